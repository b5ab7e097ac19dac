// ssu_prefill.cu -- multi-token selective state update (seq_len > 1) in one launch.
//
// Selective State Update page (TensorRT-Edge-LLM C++ API),
// mamba_ssm::invokeSelectiveStateUpdatePrefill: the decode recurrence over the tokens
// t < contextLengths[b] of a [batch, seq_len, ...] input. With the replay stash
// (replayDA, replayU, replayB, replayDT) the committed state stays read-only and the
// per-token replay inputs are written instead.
//
// The state of one (row, head) stays in registers for the whole token loop, so the pool
// is read once and (without the stash) written once; per token every state element
// costs a multiply and two FMAs, and each output row a reduction over dstate. The kernel
// is bound by FP32 issue, so the design minimises everything that is not an FMA:
//   * one CTA per (batch row, head, tile of up to 128 dim rows); a lane owns R rows x K
//     state columns (32 fp32 registers; 2 x 16 for dstate 128) in groups of 4 that
//     interleave with those of the other lanes of its row group, so a 16-byte shared load
//     of B or C serves R rows, covers consecutive addresses within the row group, and is
//     a broadcast across row groups (one wavefront per load);
//   * the update and the output partial sums use the packed two-wide FP32 instructions
//     of sm_100 (__fmul2_rn / __ffma2_rn, element-wise round-to-nearest, so each element
//     is computed exactly as by fmaf and the state matches the decode kernel bit for bit);
//   * the R partial sums of a lane are reduced across the LPR lanes sharing its rows by
//     a transposed butterfly: each step halves the values a lane holds (2 rows over 8
//     lanes take 3 shuffles);
//   * inputs are staged per chunk of TC tokens into double-buffered shared memory
//     (B and C widened to fp32, x and z, dt_eff and exp(A dt_eff)); the next chunk's raw
//     inputs are loaded into registers (as raw bits: nothing widens them before the
//     chunk ends) before the current chunk is computed, so their latency hides behind
//     TC tokens of arithmetic;
//   * per-token row sums go to shared memory, and the chunk's outputs (D skip term and
//     silu(z) gate applied) are written with coalesced stores;
//   * the replay stash is written from the staging registers (B by one CTA per group,
//     dA/dt by one CTA per head, U by every CTA for its rows);
//   * CTAs take (row, head) work in order of decreasing context length (ranked in-kernel
//     from the device lengths for batches of up to kRankMax rows, one comparison per row
//     and thread), so the longest scans start first and the tail of the launch stays
//     short; larger batches keep the natural order.
#include "ssu_common.cuh"

namespace ssu {
namespace {

constexpr int kRankMax = 32;    // batches up to this size are scheduled longest-first

// Columns of state per lane (at least N/32) and tokens per unrolled step of the scan;
// the defaults are the measured best on B200, overridable at build time for sweeps.
#ifndef SSU_PREFILL_K
#define SSU_PREFILL_K 16
#endif
#ifndef SSU_PREFILL_UNROLL
#define SSU_PREFILL_UNROLL 1
#endif
#ifndef SSU_PREFILL_PACKED
#define SSU_PREFILL_PACKED 1
#endif
constexpr int kUnroll = SSU_PREFILL_UNROLL;

template <typename S, int N> struct PGeo {
    static constexpr int KW = (N / 32) > SSU_PREFILL_K ? (N / 32) : SSU_PREFILL_K;
    static constexpr int K = KW < N ? KW : N;                // state columns per lane
    static constexpr int LPR = N / K;                        // lanes sharing a row
    static constexpr int RGW = 32 / LPR;                     // row groups per warp
    static constexpr int R = 32 / K;                         // rows per lane
    static constexpr int RPWARP = RGW * R;                   // rows per warp
    static constexpr int W = (128 / RPWARP) < 8 ? (128 / RPWARP) : 8;   // warps per CTA
    static constexpr int RTC = W * RPWARP;                   // dim rows per CTA
    static constexpr int THREADS = W * 32;
    static constexpr int TC = N > 128 ? 8 : 16;              // tokens per staged chunk
    // one staging buffer, in floats: B, C [TC][N]; x, z, row sums [TC][RTC]; dA, dt [TC]
    static constexpr int OFF_C = TC * N;
    static constexpr int OFF_X = 2 * TC * N;
    static constexpr int OFF_Z = OFF_X + TC * RTC;
    static constexpr int OFF_Y = OFF_Z + TC * RTC;
    static constexpr int OFF_DA = OFF_Y + TC * RTC;
    static constexpr int OFF_DT = OFF_DA + TC;
    static constexpr int BUF = OFF_DT + TC;
    static constexpr int SMEM = 2 * BUF * 4;
    // raw staging registers per thread: 16-byte vectors of B/C, elements of x/z
    static constexpr int VBMAX = (TC * N / 4 + THREADS - 1) / THREADS;
    static constexpr int XPT = (TC * RTC + THREADS - 1) / THREADS;
    static constexpr bool XREG = XPT <= 8;                   // else staged synchronously
    static constexpr int NVF = R >= LPR ? R / LPR : 1;       // row sums a lane ends with
    static constexpr int DUP = R >= LPR ? 1 : LPR / R;       // lanes holding the same sum
    static constexpr int XV = R % 4 == 0 ? 4 : (R % 2 == 0 ? 2 : 1);   // x floats per load
    // first column of the lane's q-th group of 4: the groups of the lanes of a row group
    // interleave, so each 16-byte shared load of B or C covers consecutive addresses
    static __device__ __forceinline__ int col(int ln, int q) { return 4 * (ln + LPR * q); }
    static_assert(K % 4 == 0 && R * K == 32 && RTC % 4 == 0 && W >= 1, "prefill geometry");
};

// Transposed butterfly over the lanes of a row group: on entry v[0..NV) are this lane's
// partial sums of NV consecutive rows; on exit v[0..) holds complete sums of the rows
// first, first+1, ... (how many: PGeo::NVF).
template <int NV, int OFF> struct Fold {
    static __device__ __forceinline__ void run(float *v, int ln, int &first)
    {
        if constexpr (OFF > 0) {
            if constexpr (NV > 1) {
                constexpr int HALF = NV / 2;
                const bool upper = (ln & OFF) != 0;
#pragma unroll
                for (int i = 0; i < HALF; ++i) {
                    const float send = upper ? v[i] : v[i + HALF];
                    const float keep = upper ? v[i + HALF] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
                }
                if (upper)
                    first += HALF;
                Fold<HALF, OFF / 2>::run(v, ln, first);
            } else {
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
                Fold<1, OFF / 2>::run(v, ln, first);
            }
        }
    }
};

__device__ __forceinline__ void widen16(const uint4 &q, int dtype, float *f)
{
    if (dtype == SSU_F32) {
        f[0] = __uint_as_float(q.x);
        f[1] = __uint_as_float(q.y);
        f[2] = __uint_as_float(q.z);
        f[3] = __uint_as_float(q.w);
    } else if (dtype == SSU_BF16) {
        Vec16<__nv_bfloat16>::unpack(q, f);
    } else {
        Vec16<__half>::unpack(q, f);
    }
}

// Length used for scheduling: padding and out-of-range rows do (almost) no work.
__device__ __forceinline__ int sched_len(const PrefillArgs &pa, int b)
{
    const int slot = pa.d.idx ? pa.d.idx[b] : b;
    if (slot < 0 || slot >= pa.d.P)
        return 0;
    const int L = pa.ctx ? pa.ctx[b] : pa.T;
    return L < 0 ? 0 : (L > pa.T ? pa.T : L);
}

template <typename S, int N>
__global__ void __launch_bounds__(PGeo<S, N>::THREADS)
ssu_prefill_kernel(const PrefillArgs pa, const int dtiles)
{
    using P = PGeo<S, N>;
    extern __shared__ __align__(16) float sm[];
    __shared__ int s_row;
    __shared__ int s_len[kRankMax];

    const DecodeArgs &a = pa.d;
    const int H = a.H, Dm = a.Dm, T = pa.T, G = a.G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---- which (row, head, dim tile): rows ranked by decreasing length
    const int per_row = H * dtiles;
    const int rank = blockIdx.x / per_row;
    const int rem = blockIdx.x % per_row;
    const int h = rem / dtiles, dtile = rem % dtiles;
    int b = rank;
    if (a.active <= kRankMax) {
        if (tid < a.active)
            s_len[tid] = sched_len(pa, tid);
        __syncthreads();
        if (tid < a.active) {
            const int mine = s_len[tid];
            int r = 0;
            for (int o = 0; o < a.active; ++o)
                r += (s_len[o] > mine) || (s_len[o] == mine && o < tid);
            if (r == rank)
                s_row = tid;
        }
        __syncthreads();
        b = s_row;
    }

    const int row0 = dtile * P::RTC;
    const bool reporter = tid == 0 && dtile == 0 && h == 0;
    const int slot = a.idx ? a.idx[b] : b;
    if (slot < 0) {                    // padding row: zero outputs at every position
        for (int i = tid; i < T * P::RTC; i += P::THREADS) {
            const int t = i / P::RTC, row = row0 + i % P::RTC;
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
    const int hpg = H / G, g = h / hpg;
    const bool write_group = stash && dtile == 0 && h % hpg == 0;
    const bool write_head = stash && dtile == 0;
    const float Ah = a.A[h];
    const float Dh = a.D ? a.D[h] : 0.f;

    // ---- this lane's rows and columns
    const int rg = lane / P::LPR, ln = lane % P::LPR;
    const int lrow = warp * P::RPWARP + rg * P::R;      // first local row of the lane
    S *base = static_cast<S *>(a.state) + (int64_t)slot * a.slot_stride + (int64_t)h * Dm * N;

    float2 st[P::R][P::K / 2];
#pragma unroll
    for (int i = 0; i < P::R; ++i) {
        const int row = row0 + lrow + i;
#pragma unroll
        for (int q = 0; q < P::K / 4; ++q) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (row < Dm)
                v = Quad<S>::load(base + (int64_t)row * N + P::col(ln, q));
            st[i][2 * q] = make_float2(v.x, v.y);
            st[i][2 * q + 1] = make_float2(v.z, v.w);
        }
    }

    // ---- staging of one chunk: raw loads into registers, then widen into a buffer
    uint4 rb[P::VBMAX], rc[P::VBMAX];
    uint32_t rx[P::XREG ? P::XPT : 1], rz[P::XREG ? P::XPT : 1];   // raw bits of x and z
    float rdt = 0.f;
    const int vb = 16 / (a.bc_dtype == SSU_F32 ? 4 : 2);   // B/C elements per 16 bytes
    const int nvec = P::TC * N / vb;

    auto load_chunk = [&](int t0) {
#pragma unroll
        for (int k = 0; k < P::VBMAX; ++k) {
            const int q = tid + k * P::THREADS;
            const int e = q * vb, t = e / N, n = e % N;
            if (q < nvec && t0 + t < L) {
                const int64_t off = (((int64_t)b * T + t0 + t) * G + g) * N + n;
                const int es = a.bc_dtype == SSU_F32 ? 4 : 2;
                rb[k] = *reinterpret_cast<const uint4 *>(static_cast<const char *>(a.B) + off * es);
                rc[k] = *reinterpret_cast<const uint4 *>(static_cast<const char *>(a.C) + off * es);
            }
        }
        if constexpr (P::XREG) {
#pragma unroll
            for (int k = 0; k < P::XPT; ++k) {
                const int e = tid + k * P::THREADS;
                const int t = e / P::RTC, row = row0 + e % P::RTC;
                rx[k] = 0u;                         // zero bits are 0.0 in every format
                rz[k] = 0u;
                if (e < P::TC * P::RTC && t0 + t < L && row < Dm) {
                    const int64_t xi = (((int64_t)b * T + t0 + t) * H + h) * Dm + row;
                    rx[k] = ld_bits(a.x, a.x_dtype, xi);
                    if (a.z)
                        rz[k] = ld_bits(a.z, a.x_dtype, xi);
                }
            }
        }
        if (tid < P::TC && t0 + tid < L)
            rdt = a.dt[((int64_t)b * T + t0 + tid) * H + h];
    };

    auto store_chunk = [&](int t0, float *buf) {
#pragma unroll
        for (int k = 0; k < P::VBMAX; ++k) {
            const int q = tid + k * P::THREADS;
            const int e = q * vb, t = e / N, n = e % N;
            if (q < nvec && t0 + t < L) {
                float fb[8], fc[8];
                widen16(rb[k], a.bc_dtype, fb);
                widen16(rc[k], a.bc_dtype, fc);
                for (int i = 0; i < vb; i += 4) {
                    const float4 b4 = make_float4(fb[i], fb[i + 1], fb[i + 2], fb[i + 3]);
                    *reinterpret_cast<float4 *>(buf + t * N + n + i) = b4;
                    *reinterpret_cast<float4 *>(buf + P::OFF_C + t * N + n + i) =
                        make_float4(fc[i], fc[i + 1], fc[i + 2], fc[i + 3]);
                    if (write_group)
                        *reinterpret_cast<float4 *>(
                            pa.st_B + (((int64_t)b * T + t0 + t) * G + g) * N + n + i) = b4;
                }
            }
        }
        for (int k = 0; k < P::XPT; ++k) {
            const int e = tid + k * P::THREADS;
            if (e >= P::TC * P::RTC)
                break;
            const int t = e / P::RTC, r = e % P::RTC, row = row0 + r;
            float xv = 0.f, zv = 0.f;
            const bool in = t0 + t < L && row < Dm;
            const int64_t xi = (((int64_t)b * T + t0 + t) * H + h) * Dm + row;
            if constexpr (P::XREG) {
                xv = bits_f32(rx[k], a.x_dtype);
                zv = bits_f32(rz[k], a.x_dtype);
            } else if (in) {
                xv = ld_f32(a.x, a.x_dtype, xi);
                if (a.z)
                    zv = ld_f32(a.z, a.x_dtype, xi);
            }
            buf[P::OFF_X + t * P::RTC + r] = xv;
            buf[P::OFF_Z + t * P::RTC + r] = zv;
            if (stash && in)
                pa.st_U[xi] = xv;
        }
        if (tid < P::TC && t0 + tid < L) {
            const int64_t bth = ((int64_t)b * T + t0 + tid) * H + h;
            const float dte = effective_dt(rdt, a.dt_bias, h, a.softplus);
            const float dA = expf(Ah * dte);
            buf[P::OFF_DT + tid] = dte;
            buf[P::OFF_DA + tid] = dA;
            if (write_head) {
                pa.st_dA[bth] = dA;
                pa.st_dt[bth] = dte;
            }
        }
    };

    load_chunk(0);
    store_chunk(0, sm);
    __syncthreads();

    for (int c = 0, t0 = 0; t0 < L; ++c, t0 += P::TC) {
        float *cur = sm + (c & 1) * P::BUF;
        float *nxt = sm + ((c & 1) ^ 1) * P::BUF;
        const int nt = min(P::TC, L - t0);
        const bool more = t0 + P::TC < L;
        if (more)
            load_chunk(t0 + P::TC);            // in flight during this chunk's arithmetic

        // ---- the recurrence, token by token, state in registers
        auto token = [&](const int t) {
            const float dA = cur[P::OFF_DA + t];
            const float dte = cur[P::OFF_DT + t];
            const float2 dA2 = make_float2(dA, dA);
            float2 B2[P::K / 2], C2[P::K / 2];
#pragma unroll
            for (int q = 0; q < P::K / 4; ++q) {
                const float4 b4 = *reinterpret_cast<const float4 *>(cur + t * N + P::col(ln, q));
                const float4 c4 =
                    *reinterpret_cast<const float4 *>(cur + P::OFF_C + t * N + P::col(ln, q));
                B2[2 * q] = make_float2(b4.x, b4.y);
                B2[2 * q + 1] = make_float2(b4.z, b4.w);
                C2[2 * q] = make_float2(c4.x, c4.y);
                C2[2 * q + 1] = make_float2(c4.z, c4.w);
            }
            float xv[P::R];
            const float *xt = cur + P::OFF_X + t * P::RTC + lrow;
#pragma unroll
            for (int q = 0; q < P::R; q += P::XV) {
                if constexpr (P::XV == 4) {
                    const float4 x4 = *reinterpret_cast<const float4 *>(xt + q);
                    xv[q] = x4.x;
                    xv[q + 1] = x4.y;
                    xv[q + 2] = x4.z;
                    xv[q + 3] = x4.w;
                } else if constexpr (P::XV == 2) {
                    const float2 x2 = *reinterpret_cast<const float2 *>(xt + q);
                    xv[q] = x2.x;
                    xv[q + 1] = x2.y;
                } else {
                    xv[q] = xt[q];
                }
            }
            float part[P::R];
#pragma unroll
            for (int i = 0; i < P::R; ++i) {
                const float dtx = dte * xv[i];
                const float2 d2 = make_float2(dtx, dtx);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < P::K / 2; ++k) {
#if SSU_PREFILL_PACKED
                    st[i][k] = __ffma2_rn(st[i][k], dA2, __fmul2_rn(B2[k], d2));
                    acc = __ffma2_rn(st[i][k], C2[k], acc);
#else
                    st[i][k].x = fmaf(st[i][k].x, dA, B2[k].x * dtx);
                    st[i][k].y = fmaf(st[i][k].y, dA, B2[k].y * dtx);
                    acc.x = fmaf(st[i][k].x, C2[k].x, acc.x);
                    acc.y = fmaf(st[i][k].y, C2[k].y, acc.y);
#endif
                }
                part[i] = acc.x + acc.y;
            }
            int first = 0;
            Fold<P::R, P::LPR / 2>::run(part, ln, first);
            if (ln % P::DUP == 0) {
#pragma unroll
                for (int i = 0; i < P::NVF; ++i)
                    cur[P::OFF_Y + t * P::RTC + lrow + first + i] = part[i];
            }
        };
        int t = 0;
        for (; t + kUnroll <= nt; t += kUnroll) {
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                token(t + u);
        }
        for (; t < nt; ++t)
            token(t);
        __syncthreads();                         // row sums of this chunk complete

        // ---- outputs of the chunk: skip term and gate, coalesced along dim
        for (int i = tid; i < nt * P::RTC; i += P::THREADS) {
            const int t = i / P::RTC, r = i % P::RTC, row = row0 + r;
            if (row < Dm) {
                float y = cur[P::OFF_Y + t * P::RTC + r] + Dh * cur[P::OFF_X + t * P::RTC + r];
                if (a.z)
                    y *= silu_f(cur[P::OFF_Z + t * P::RTC + r]);
                st_f32(a.out, a.x_dtype, (((int64_t)b * T + t0 + t) * H + h) * Dm + row, y);
            }
        }
        if (more)
            store_chunk(t0 + P::TC, nxt);
        __syncthreads();                         // next chunk staged; this one consumed
    }

    // ---- final state, once (the stash mode leaves the committed state read-only)
    if (!stash) {
#pragma unroll
        for (int i = 0; i < P::R; ++i) {
            const int row = row0 + lrow + i;
            if (row < Dm) {
#pragma unroll
                for (int q = 0; q < P::K / 4; ++q)
                    Quad<S>::store(base + (int64_t)row * N + P::col(ln, q),
                                   make_float4(st[i][2 * q].x, st[i][2 * q].y,
                                               st[i][2 * q + 1].x, st[i][2 * q + 1].y));
            }
        }
    }
}

template <typename S, int N>
int launch_n(const PrefillArgs &a, cudaStream_t s)
{
    using P = PGeo<S, N>;
    const int64_t dtiles = (a.d.Dm + P::RTC - 1) / P::RTC;
    const int64_t grid = (int64_t)a.d.active * a.d.H * dtiles;
    if (grid == 0 || a.T == 0)
        return SSU_OK;
    if (grid > 0x7fffffffLL)
        return SSU_ERR_SHAPE;
    static bool configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        dev = 0;
    if (!configured[dev]) {
        cudaFuncSetAttribute(ssu_prefill_kernel<S, N>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM);
        configured[dev] = true;
    }
    ssu_prefill_kernel<S, N><<<(unsigned)grid, P::THREADS, P::SMEM, s>>>(a, (int)dtiles);
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
