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
// costs a multiply and two FMAs. The kernel is bound by FP32 issue, so the design spends
// as few instructions as possible on anything else:
//   * a lane owns whole state rows (all N columns of R rows, 128 fp32 registers at
//     dstate 128; above 128 columns two lanes share a row). The dstate reduction of an
//     output row then completes inside the lane -- no shuffles -- and every lane of a
//     warp reads the same B and C values, so each 16-byte shared load is a broadcast
//     (one wavefront);
//   * the update and the output sums use the packed two-wide FP32 instructions of sm_100
//     (__fmul2_rn / __ffma2_rn, element-wise round-to-nearest, so every element is
//     computed exactly as fmaf(s, dA, B * (dt * x)) and the state matches the decode
//     kernel bit for bit), with four partial sums per row to shorten dependency chains;
//   * inputs arrive per chunk of kTC tokens: B, C, x and z are fetched by the bulk-copy
//     engine (cp.async.bulk, completion on an mbarrier, bounded waits) into a
//     double-buffered raw stage one chunk ahead; B and C are widened to fp32 once per
//     chunk; x and z are widened where they are used; shapes whose rows are not 16-byte
//     aligned take a plain-load path instead;
//   * outputs (D skip term and silu(z) gate applied) and the U stash are written by the
//     lane that owns the row, 32 consecutive rows per warp store;
//   * CTAs of two warps with a register budget that keeps several CTAs per SM resident,
//     so each scheduler has more than one warp of FMAs to interleave;
//   * CTAs take (row, head) work in order of decreasing context length (ranked in-kernel
//     from the device lengths for batches of up to kRankMax rows), so the longest scans
//     start first.
#include "ssu_async.cuh"
#include "ssu_common.cuh"

namespace ssu {
namespace {

// Tokens per staged chunk and the register budget (CTAs of kWarpsPerCta warps that must
// fit kMinCtas per SM); the defaults are the measured best on B200, overridable at build
// time for tuning sweeps.
#ifndef SSU_PREFILL_TC
#define SSU_PREFILL_TC 16
#endif
#ifndef SSU_PREFILL_MIN_CTAS
#define SSU_PREFILL_MIN_CTAS 4
#endif
#ifndef SSU_PREFILL_NA
#define SSU_PREFILL_NA 4
#endif
#ifndef SSU_PREFILL_UNROLL_T
#define SSU_PREFILL_UNROLL_T 1
#endif
#define SSU_STRINGIFY(x) #x
#define SSU_PRAGMA_UNROLL(n) _Pragma(SSU_STRINGIFY(unroll n))
constexpr int kTC = SSU_PREFILL_TC;
constexpr int kWarpsPerCta = 2;
constexpr int kMinCtas = SSU_PREFILL_MIN_CTAS;

template <int N> struct PGeo {
    static constexpr int LPR = N > 128 ? N / 128 : 1;        // lanes sharing a row
    static constexpr int K = N / LPR;                        // state columns per lane
    static constexpr int R = N >= 128 ? 1 : ((128 / N) < 4 ? (128 / N) : 4);   // rows/lane
    static constexpr int RSTEP = 32 / LPR;                   // row stride inside a warp
    static constexpr int RW = RSTEP * R;                     // rows per warp
    static constexpr int NA = SSU_PREFILL_NA < K / 4 ? SSU_PREFILL_NA : K / 4;  // partial sums
    static_assert(K % 4 == 0 && (K / 4) % NA == 0, "prefill geometry");
};

// Shared-memory layout of one CTA, all offsets 16-byte aligned: two raw stages (B, C, x,
// z in their storage types), B and C widened to fp32, dA and dt_eff per token, barriers.
struct PLayout {
    int raw_b, raw_c, raw_x, raw_z, raw_bytes;
    int f_b, f_c, f_da, f_dt, bars, total;
    __host__ __device__ static int up16(int v) { return (v + 15) & ~15; }
    __host__ __device__ PLayout(int N, int rtc, int es_bc, int es_x)
    {
        raw_b = 0;
        raw_c = up16(kTC * N * es_bc);
        raw_x = raw_c + up16(kTC * N * es_bc);
        raw_z = raw_x + up16(kTC * rtc * es_x);
        raw_bytes = raw_z + up16(kTC * rtc * es_x);
        f_b = 2 * raw_bytes;
        f_c = f_b + kTC * N * 4;
        f_da = f_c + kTC * N * 4;
        f_dt = f_da + kTC * 4;
        bars = up16(f_dt + kTC * 4);
        total = bars + 16;
    }
};

template <typename S, int N>
__global__ void __launch_bounds__(kWarpsPerCta * 32, kMinCtas)
ssu_prefill_kernel(const PrefillArgs pa, const int dtiles, const int rtc, const int bulk)
{
    using P = PGeo<N>;
    extern __shared__ __align__(16) uint8_t sm[];
    __shared__ int s_row;
    __shared__ int s_len[kRankMax];

    const DecodeArgs &a = pa.d;
    const int H = a.H, Dm = a.Dm, T = pa.T, G = a.G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthreads = blockDim.x;
    const int es_bc = a.bc_dtype == SSU_F32 ? 4 : 2;
    const int es_x = a.x_dtype == SSU_F32 ? 4 : 2;
    const PLayout lay(N, rtc, es_bc, es_x);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + lay.bars);
    float *fB = reinterpret_cast<float *>(sm + lay.f_b);
    float *fC = reinterpret_cast<float *>(sm + lay.f_c);
    float *sdA = reinterpret_cast<float *>(sm + lay.f_da);
    float *sdt = reinterpret_cast<float *>(sm + lay.f_dt);

    // ---- which (row, head, dim tile): rows ranked by decreasing length
    const int per_row = H * dtiles;
    const int rank = blockIdx.x / per_row;
    const int rem = blockIdx.x % per_row;
    const int h = rem / dtiles, dtile = rem % dtiles;
    const int b = prefill_ranked_row(pa, rank, s_len, &s_row);

    const int row0 = dtile * rtc;
    const int rows_c = min(rtc, Dm - row0);
    const bool reporter = tid == 0 && dtile == 0 && h == 0;
    const int slot = a.idx ? a.idx[b] : b;
    if (slot < 0) {                    // padding row: zero outputs at every position
        for (int i = tid; i < T * rows_c; i += nthreads) {
            const int t = i / rows_c, row = row0 + i % rows_c;
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
    const char *Bg = static_cast<const char *>(a.B);
    const char *Cg = static_cast<const char *>(a.C);
    const char *Xg = static_cast<const char *>(a.x);
    const char *Zg = static_cast<const char *>(a.z);

    // ---- fetch chunk c (tokens c*kTC ..) into raw stage c & 1
    auto fetch = [&](int c) {
        uint8_t *raw = sm + (c & 1) * lay.raw_bytes;
        const int t0 = c * kTC, nt = min(kTC, L - t0);
        const int64_t bt0 = (int64_t)b * T + t0;
        if (bulk) {                    // one thread drives the copy engine
            if (tid == 0) {
                uint64_t *bar = &full[c & 1];
                const uint32_t nb = (uint32_t)(N * es_bc), nx = (uint32_t)(rows_c * es_x);
                mbar_arrive_expect_tx(bar, 2u * nt * nb + (a.z ? 2u : 1u) * nt * nx +
                                               fault_tx(kFaultPrefill, -1, c));
                if (G == 1) {
                    bulk_load(raw + lay.raw_b, Bg + bt0 * nb, nt * nb, bar);
                    bulk_load(raw + lay.raw_c, Cg + bt0 * nb, nt * nb, bar);
                } else {
                    for (int t = 0; t < nt; ++t) {
                        const int64_t off = ((bt0 + t) * G + g) * nb;
                        bulk_load(raw + lay.raw_b + t * nb, Bg + off, nb, bar);
                        bulk_load(raw + lay.raw_c + t * nb, Cg + off, nb, bar);
                    }
                }
                for (int t = 0; t < nt; ++t) {
                    const int64_t off = (((bt0 + t) * H + h) * Dm + row0) * es_x;
                    bulk_load(raw + lay.raw_x + t * rtc * es_x, Xg + off, nx, bar);
                    if (a.z)
                        bulk_load(raw + lay.raw_z + t * rtc * es_x, Zg + off, nx, bar);
                }
            }
        } else {                       // rows not 16-byte aligned: plain loads, synchronous
            for (int i = tid; i < nt * N; i += nthreads) {
                const int t = i / N, n = i % N;
                const int64_t off = ((bt0 + t) * G + g) * N + n;
                memcpy(raw + lay.raw_b + (t * N + n) * es_bc, Bg + off * es_bc, es_bc);
                memcpy(raw + lay.raw_c + (t * N + n) * es_bc, Cg + off * es_bc, es_bc);
            }
            for (int i = tid; i < nt * rows_c; i += nthreads) {
                const int t = i / rows_c, r = i % rows_c;
                const int64_t off = ((bt0 + t) * H + h) * Dm + row0 + r;
                memcpy(raw + lay.raw_x + (t * rtc + r) * es_x, Xg + off * es_x, es_x);
                if (a.z)
                    memcpy(raw + lay.raw_z + (t * rtc + r) * es_x, Zg + off * es_x, es_x);
            }
        }
    };

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        fence_mbar_init();
    }
    __syncthreads();

    // ---- this lane's rows and columns: rows rbase + i*RSTEP, float4 groups q*LPR + ln
    const int ln = lane % P::LPR;
    const int rbase = warp * P::RW + lane / P::LPR;
    S *base = static_cast<S *>(a.state) + (int64_t)slot * a.slot_stride + (int64_t)h * Dm * N;
    float2 st[P::R][P::K / 2];
#pragma unroll
    for (int i = 0; i < P::R; ++i) {
        const int r = rbase + i * P::RSTEP;
        const bool in = r < rows_c;
#pragma unroll
        for (int q = 0; q < P::K / 4; ++q) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (in)
                v = Quad<S>::load(base + (int64_t)(row0 + r) * N + 4 * (q * P::LPR + ln));
            st[i][2 * q] = make_float2(v.x, v.y);
            st[i][2 * q + 1] = make_float2(v.z, v.w);
        }
    }

    const int nchunks = (L + kTC - 1) / kTC;
    fetch(0);
    if (nchunks > 1)
        fetch(1);
    float rdt = 0.f;                                     // dt of the coming chunk (tid < kTC)
    if (tid < kTC && tid < L)
        rdt = a.dt[((int64_t)b * T + tid) * H + h];
    const int ve = 16 / es_bc;                           // B/C elements per 16 bytes

    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * kTC, nt = min(kTC, L - t0);
        const uint8_t *raw = sm + (c & 1) * lay.raw_bytes;
        if (bulk) {
            if (!__syncthreads_and(mbar_wait(&full[c & 1], (uint32_t)(c >> 1) & 1u))) {
                // Never expected: report, wait (bounded) for both chunks in flight so
                // that their copies land before the CTA ends, stop.
                if (tid == 0) {
                    if (a.err)
                        atomicOr(a.err, SSU_FLAG_TIMEOUT);
                    for (int cc = c; cc < min(c + 2, nchunks); ++cc)
                        mbar_wait(&full[cc & 1], (uint32_t)(cc >> 1) & 1u);
                }
                return;
            }
        } else {
            __syncthreads();
        }
        // ---- widen B and C (16 bytes at a time), finish dt and dA, write the token stash
        for (int i = tid * ve; i < nt * N; i += nthreads * ve) {
            float fb[8], fc[8];
            const uint4 qb = *reinterpret_cast<const uint4 *>(raw + lay.raw_b + i * es_bc);
            const uint4 qc = *reinterpret_cast<const uint4 *>(raw + lay.raw_c + i * es_bc);
            if (a.bc_dtype == SSU_F32) {
                Vec16<float>::unpack(qb, fb);
                Vec16<float>::unpack(qc, fc);
            } else if (a.bc_dtype == SSU_BF16) {
                Vec16<__nv_bfloat16>::unpack(qb, fb);
                Vec16<__nv_bfloat16>::unpack(qc, fc);
            } else {
                Vec16<__half>::unpack(qb, fb);
                Vec16<__half>::unpack(qc, fc);
            }
            for (int e = 0; e < ve; e += 4) {
                const float4 b4 = make_float4(fb[e], fb[e + 1], fb[e + 2], fb[e + 3]);
                *reinterpret_cast<float4 *>(fB + i + e) = b4;
                *reinterpret_cast<float4 *>(fC + i + e) =
                    make_float4(fc[e], fc[e + 1], fc[e + 2], fc[e + 3]);
                if (write_group)
                    *reinterpret_cast<float4 *>(
                        pa.st_B + (((int64_t)b * T + t0 + (i + e) / N) * G + g) * N +
                        (i + e) % N) = b4;
            }
        }
        if (tid < nt) {
            const int64_t bth = ((int64_t)b * T + t0 + tid) * H + h;
            const float dte = effective_dt(rdt, a.dt_bias, h, a.softplus);
            const float dA = expf(Ah * dte);
            sdt[tid] = dte;
            sdA[tid] = dA;
            if (write_head) {
                pa.st_dA[bth] = dA;
                pa.st_dt[bth] = dte;
            }
            if (t0 + kTC + tid < L)                      // prefetch the next chunk's dt
                rdt = a.dt[((int64_t)b * T + t0 + kTC + tid) * H + h];
        }
        __syncthreads();

        // ---- the recurrence, token by token, state in registers
        SSU_PRAGMA_UNROLL(SSU_PREFILL_UNROLL_T)
        for (int t = 0; t < nt; ++t) {
            const float dA = sdA[t];
            const float dte = sdt[t];
            const float2 dA2 = make_float2(dA, dA);
            float xv[P::R];
            float2 d2[P::R];
            float2 acc[P::R][P::NA];
#pragma unroll
            for (int i = 0; i < P::R; ++i) {
                const int r = rbase + i * P::RSTEP;
                xv[i] = r < rows_c ? ld_f32(raw + lay.raw_x, a.x_dtype, t * rtc + r) : 0.f;
                const float dtx = dte * xv[i];
                d2[i] = make_float2(dtx, dtx);
#pragma unroll
                for (int j = 0; j < P::NA; ++j)
                    acc[i][j] = make_float2(0.f, 0.f);
            }
            const float *Bt = fB + t * N;
            const float *Ct = fC + t * N;
#pragma unroll
            for (int q = 0; q < P::K / 4; ++q) {
                const float4 b4 = *reinterpret_cast<const float4 *>(Bt + 4 * (q * P::LPR + ln));
                const float4 c4 = *reinterpret_cast<const float4 *>(Ct + 4 * (q * P::LPR + ln));
                const float2 b01 = make_float2(b4.x, b4.y), b23 = make_float2(b4.z, b4.w);
                const float2 c01 = make_float2(c4.x, c4.y), c23 = make_float2(c4.z, c4.w);
#pragma unroll
                for (int i = 0; i < P::R; ++i) {
                    st[i][2 * q] = __ffma2_rn(st[i][2 * q], dA2, __fmul2_rn(b01, d2[i]));
                    st[i][2 * q + 1] = __ffma2_rn(st[i][2 * q + 1], dA2, __fmul2_rn(b23, d2[i]));
                    acc[i][q % P::NA] = __ffma2_rn(st[i][2 * q], c01, acc[i][q % P::NA]);
                    acc[i][q % P::NA] = __ffma2_rn(st[i][2 * q + 1], c23, acc[i][q % P::NA]);
                }
            }
#pragma unroll
            for (int i = 0; i < P::R; ++i) {
                float y = 0.f;
#pragma unroll
                for (int j = 0; j < P::NA; ++j)
                    y += acc[i][j].x + acc[i][j].y;
                if constexpr (P::LPR > 1)
                    y += __shfl_xor_sync(0xffffffffu, y, 1);
                const int r = rbase + i * P::RSTEP;
                if (ln == 0 && r < rows_c) {
                    const int64_t xi = (((int64_t)b * T + t0 + t) * H + h) * Dm + row0 + r;
                    y += Dh * xv[i];
                    if (a.z) {
                        // silu(z) = z * sigmoid(z), with the fast exponential and division
                        // (relative error ~1e-7, far inside the output tolerance)
                        const float zv = ld_f32(raw + lay.raw_z, a.x_dtype, t * rtc + r);
                        y *= __fdividef(zv, 1.f + __expf(-zv));
                    }
                    st_f32(a.out, a.x_dtype, xi, y);
                    if (stash)
                        pa.st_U[xi] = xv[i];
                }
            }
        }
        __syncthreads();                                 // raw stage c & 1 and fB/fC free
        if (c + 2 < nchunks)
            fetch(c + 2);
    }

    // ---- final state, once (the stash mode leaves the committed state read-only)
    if (!stash) {
#pragma unroll
        for (int i = 0; i < P::R; ++i) {
            const int r = rbase + i * P::RSTEP;
            if (r < rows_c) {
#pragma unroll
                for (int q = 0; q < P::K / 4; ++q)
                    Quad<S>::store(base + (int64_t)(row0 + r) * N + 4 * (q * P::LPR + ln),
                                   make_float4(st[i][2 * q].x, st[i][2 * q].y,
                                               st[i][2 * q + 1].x, st[i][2 * q + 1].y));
            }
        }
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Shared memory of the largest prefill layout at dstate N (fp32 B/C, x and z).
template <int N>
int smem_limit()
{
    return PLayout(N, kWarpsPerCta * PGeo<N>::RW, 4, 4).total;
}

template <typename S, int N>
int launch_n(const PrefillArgs &a, cudaStream_t s)
{
    using P = PGeo<N>;
    const int Dm = a.d.Dm;
    const int warps = kWarpsPerCta;
    const int rtc = warps * P::RW;
    const int64_t dtiles = (Dm + rtc - 1) / rtc;
    const int64_t grid = (int64_t)a.d.active * a.d.H * dtiles;
    if (grid == 0 || a.T == 0)
        return SSU_OK;
    if (grid > 0x7fffffffLL)
        return SSU_ERR_SHAPE;
    const int es_bc = a.d.bc_dtype == SSU_F32 ? 4 : 2;
    const int es_x = a.d.x_dtype == SSU_F32 ? 4 : 2;
    // Bulk copies need 16-byte aligned rows: B/C rows always are (N >= 8 elements of at
    // least 2 bytes, 16-byte aligned base checked by the caller); x/z rows are when Dm
    // and the dim tile are multiples of 16 bytes.
    const int bulk = aligned16(a.d.x) && (!a.d.z || aligned16(a.d.z)) &&
                     (Dm * es_x) % 16 == 0 && (rtc * es_x) % 16 == 0;
    const PLayout lay(N, rtc, es_bc, es_x);
    // the limit is raised once to the largest layout any dtype combination needs
    const KernelFacts *f = kernel_facts<ssu_prefill_kernel<S, N>>(warps * 32, smem_limit<N>());
    if (!f || f->status != SSU_OK || lay.total > smem_limit<N>())
        return SSU_ERR_CUDA;
    return launch_kernel(ssu_prefill_kernel<S, N>, (unsigned)grid, warps * 32, lay.total, s, a,
                         (int)dtiles, rtc, bulk);
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

#ifdef SSU_WAIT_TEST
SSU_WAIT_FAULT_SETTER(wait_fault_set_prefill)
#endif

int launch_prefill(const PrefillArgs &a, int state_dtype, cudaStream_t s)
{
    const int tc = launch_prefill_tc(a, state_dtype, s);   // the chunked tensor-core form
    if (tc >= 0)
        return tc;
    switch (state_dtype) {
    case SSU_F32: return launch_s<float>(a, s);
    case SSU_F16: return launch_s<__half>(a, s);
    case SSU_BF16: return launch_s<__nv_bfloat16>(a, s);
    default: return SSU_ERR_DTYPE;
    }
}

}  // namespace ssu
