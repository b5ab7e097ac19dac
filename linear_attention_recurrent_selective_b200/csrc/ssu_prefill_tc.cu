// ssu_prefill_tc.cu -- the multi-token prefill on the tcgen05 tensor cores (chunked form).
//
// Selective State Update page (TensorRT-Edge-LLM C++ API),
// mamba_ssm::invokeSelectiveStateUpdatePrefill: the decode recurrence
//     s_t = a_t s_{t-1} + dt_t x_t B_t^T,   y_t = s_t C_t + D x_t  (times silu(z_t)),
//     a_t = exp(A dt_t),
// over the tokens t < contextLengths[b] of one launch, with the optional replay stash. The
// contract is the one of ssu_prefill.cu; this file evaluates the same recurrence in another
// order. Over a chunk of up to L = 128 tokens, with Lambda_t = sum over l <= t of A dt_l
// (counted from the chunk's start, in double) and w(t, m) = exp(Lambda_t - Lambda_m), the
// product of the decays of tokens m+1 .. t, the state s at the chunk's start unrolls to
//     y_t   = e^{Lambda_t} (C_t . s) + sum_{m <= t} w(t, m) dt_m (C_t . B_m) x_m + D x_t
//     s_end = e^{Lambda_last} s + sum_m w(last, m) dt_m x_m B_m^T
// whose dense parts are four matrix products per (row, head, 64-row dim tile) and chunk,
// each a chain of tcgen05.mma (kind::f16, bf16 operands from shared memory in the
// K-major 128-byte-swizzled layout, fp32 accumulators in tensor memory):
//     D1[t][d] = sum_n C[t][n] s[d][n]              A = C, B = s in three bf16 pieces
//     D2[t][m] = sum_n C[t][n] B[m][n]              A = C, B = B
//     D3[t][d] = sum_m G[t][m] X[m][d]              A = G in three bf16 pieces, B = X^T
//         with G[t][m] = D2[t][m] w(t, m) dt_m for m <= t, else 0
//     D4[n][d] = sum_m B[m][n] w(last, m) dt_m X[m][d]   A = B^T, B = (w dt X)^T in pieces
// after which y = e^{Lambda_t} D1 + D3 + D x (gated) and s_end = e^{Lambda_last} s + D4^T.
// Every fp32 operand (the state, G, w dt X) is split into three bf16 pieces that sum to it
// exactly (p1 = v with its low 16 bits cleared, p2 the same of v - p1, p3 = v - p1 - p2:
// each difference exact in fp32, p3 within the 8 significant bits of a bf16); bf16 inputs
// enter exactly; products of two bf16 values are exact in the fp32 accumulator. Where the
// pieces are the B operand (D1, D4) they are stacked as one operand of 192 rows, so one
// chain of N = 192 gives the three partial products side by side; G's pieces, the A
// operand of D3, take a chain each. The results therefore carry fp32 accuracy: the same
// values as the sequential form up to the order of the fp32 sums. (Two pieces, 2^-17, were
// measured not to be enough even for the bf16 outputs: the error is relative to the terms
// summed, and where terms of order 10 cancel to an output near zero it exceeds the 1e-5
// absolute part of the tolerance.)
//
// Work: one CTA of 8 warps per (row, head, dim tile), rows ranked longest first; the
// state lives in registers (thread (n, half) holds s[d][n] for 32 dim rows d) and in
// shared memory as the three pieces of the next D1. Per chunk: the chunk's C, B and x rows
// arrive by cp.async (issued while the previous chunk's epilogue runs); one thread issues
// D1 and D2 while the others transpose B and x into B^T and X^T; G and (w dt X)^T are
// formed over the buffers the first products no longer need; one thread issues D3 and D4;
// then every thread finishes its token's outputs and its state column. Shared memory is
// reused across the phases (C and B, then G; the state pieces, then (w dt X)^T), 211 KB
// in all, one CTA per SM holding the whole tensor memory.
//
// Applies to bf16 x (and z), bf16 B and C, dstate 128 and dim a multiple of 8 with
// 16-byte aligned rows; every other case runs the CUDA-core form of ssu_prefill.cu.
#include "ssu_async.cuh"
#include "ssu_common.cuh"
#include "ssu_tc.cuh"

namespace ssu {
namespace {

constexpr int kL = 128;                 // tokens per chunk: M of every product
constexpr int kDT = 64;                 // dim rows per CTA: N of D1, D3, D4
constexpr int kNS = 128;                // dstate
constexpr int kThr = 256;               // 8 warps; warp w reads TMEM lanes 32 (w % 4) ..
constexpr uint32_t kCols = 512;         // tensor-memory columns, the whole SM's
// Accumulator columns. D1 and D4 take the three pieces of their B operand stacked as one
// operand of 192 rows (64 per piece), so each is one MMA chain of N = 192 whose three
// 64-column blocks are summed in the epilogue; D4 reuses D2's columns, which phase 2 has
// read before phase 3 issues it.
constexpr uint32_t kD1 = 0, kD3 = 192, kD2 = 256, kD4 = 256;

// bf16 pieces per operand (G, the state's copy in D1, (w dt X)^T)
constexpr int kPG = 3, kPS = 3, kPW = 3;

// Shared memory, byte offsets from a 1024-byte aligned base. A K-block (64 columns) of a
// 128-row bf16 operand is kBlkM bytes, of a 64-row one kBlkN.
constexpr int kBlkM = kL * 128;
constexpr int kBlkN = kDT * 128;
constexpr int kOffC = 0;                          // C chunk [t][n]            (phase 1)
constexpr int kOffB = kOffC + 2 * kBlkM;          // B chunk [m][n]            (phase 1)
constexpr int kOffG = 0;                          // G pieces [t][m]           (phase 2)
constexpr int kPieceG = 2 * kBlkM;
constexpr int kOffS = kOffG + kPG * kPieceG;      // state pieces [d][n]       (phase 1)
constexpr int kOffW = kOffS;                      // (w dt X)^T pieces [d][m]  (phase 2)
constexpr int kPieceN = 2 * kBlkN;
constexpr int kOffBT = kOffS + kPW * kPieceN;     // B^T [n][m]
constexpr int kOffXT = kOffBT + 2 * kBlkM;        // X^T [d][m]
constexpr int kOffX = kOffXT + kPieceN;           // x rows [t][d], 128 B a row (epilogue;
                                                   // chunks swizzled by t % 8)
constexpr int kOffXL = kOffG + 2 * kPieceG;       // where the next chunk's x rows land: in
                                                  // the third G piece, free from the last
                                                  // products' completion to phase 2
constexpr int kOffLam = kOffX + kL * kDT * 2;     // Lambda_t (log2 units) as a float pair
constexpr int kOffDt = kOffLam + kL * 8;          // dt_eff of each token
constexpr int kOffPt = kOffDt + kL * 4;           // e^{Lambda_t}
constexpr int kOffWl = kOffPt + kL * 4;           // w(last, m) dt_m
constexpr int kOffTot = kOffWl + kL * 4;          // per-warp Lambda totals (4 doubles)
static_assert(kPG * kPieceG >= kOffB + 2 * kBlkM && kPS <= kPW, "G over C and B");
constexpr int kOffBar = kOffTot + 32;             // two mbarriers: D1 and D2, D3 and D4
constexpr int kOffTptr = kOffBar + 16;
constexpr int kSmem = kOffTptr + 16 + 1024;       // + slack for aligning the base
constexpr double kLog2e = 1.4426950408889634;
static_assert(kOffS % 1024 == 0 && kOffBT % 1024 == 0 && kOffXT % 1024 == 0,
              "operands start on 1024-byte boundaries");
static_assert(kSmem <= 227 * 1024, "shared memory of the chunked prefill");

__device__ __forceinline__ void zero16(uint8_t *p)
{
    *reinterpret_cast<uint4 *>(p) = make_uint4(0u, 0u, 0u, 0u);
}

// 8 x 8 transpose of 16-bit values: in[i] is row i (8 values), out[j] is column j.
__device__ __forceinline__ void transpose8(const uint4 (&in)[8], uint4 (&out)[8])
{
    uint32_t a[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        a[i][0] = in[i].x;
        a[i][1] = in[i].y;
        a[i][2] = in[i].z;
        a[i][3] = in[i].w;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t o[4];
#pragma unroll
        for (int w = 0; w < 4; ++w)
            o[w] = __byte_perm(a[2 * w][j >> 1], a[2 * w + 1][j >> 1],
                               (j & 1) ? 0x7632 : 0x5410);
        out[j] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// NP bf16 pieces of eight fp32 values, packed 16 bytes each. Each piece is the rest so
// far with its low 16 bits cleared (bf16 truncation), and the rest after it is exact (the
// cleared bits); three pieces hold an fp32 value exactly.
template <int NP>
__device__ __forceinline__ void split8(const float (&v)[8], uint4 (&p)[NP])
{
    float r[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        r[e] = v[e];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t u0 = __float_as_uint(r[2 * q]), u1 = __float_as_uint(r[2 * q + 1]);
            w[q] = __byte_perm(u0, u1, 0x7632);      // the two high halves
            if (k + 1 < NP) {
                r[2 * q] -= __uint_as_float(u0 & 0xFFFF0000u);
                r[2 * q + 1] -= __uint_as_float(u1 & 0xFFFF0000u);
            }
        }
        p[k] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// 2^v by the special-function unit (ex2.approx.ftz: about 2^-22 relative error, results
// below 2^-126 flushed to zero, which is what a decay that small contributes anyway).
__device__ __forceinline__ float pow2(float v)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

// The ssu_dtype code of a state storage type.
template <typename S> struct StateCode { static constexpr int v = SSU_F32; };
template <> struct StateCode<__half> { static constexpr int v = SSU_F16; };
template <> struct StateCode<__nv_bfloat16> { static constexpr int v = SSU_BF16; };

// NP bf16 pieces of one fp32 value (truncation, as split8).
template <int NP>
__device__ __forceinline__ void split1(float v, __nv_bfloat16 (&p)[NP])
{
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const uint32_t u = __float_as_uint(v);
        p[k] = __ushort_as_bfloat16(static_cast<unsigned short>(u >> 16));
        v -= __uint_as_float(u & 0xFFFF0000u);
    }
}

template <typename S>
__global__ void __launch_bounds__(kThr, 1)
ssu_prefill_tc_kernel(const __grid_constant__ PrefillArgs pa, const int dtiles)
{
    extern __shared__ __align__(16) uint8_t sm_dyn[];
    uint8_t *sm = sm_dyn + ((1024 - (smem_u32(sm_dyn) & 1023)) & 1023);
    __shared__ int s_row;
    __shared__ int s_len[kRankMax];

    const DecodeArgs &a = pa.d;
    const int H = a.H, Dm = a.Dm, T = pa.T, G = a.G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, half = warp >> 2;
    const int r = 32 * quarter + lane;    // this thread's TMEM lane: token t, or state column n

    // ---- which (row, head, dim tile)
    const int per_row = H * dtiles;
    const int rank = blockIdx.x / per_row;
    const int h = (blockIdx.x % per_row) / dtiles, dtile = blockIdx.x % dtiles;
    const int b = prefill_ranked_row(pa, rank, s_len, &s_row);
    const int row0 = dtile * kDT, rows = min(kDT, Dm - row0);
    const bool reporter = tid == 0 && dtile == 0 && h == 0;
    const int slot = a.idx ? a.idx[b] : b;
    if (slot < 0) {                          // padding row: zero outputs at every position
        for (int i = tid; i < T * rows; i += kThr) {
            const int t = i / rows, d = row0 + i % rows;
            st_f32(a.out, a.x_dtype, (((int64_t)b * T + t) * H + h) * Dm + d, 0.f);
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
    const __nv_bfloat16 *Cg = static_cast<const __nv_bfloat16 *>(a.C);
    const __nv_bfloat16 *Bg = static_cast<const __nv_bfloat16 *>(a.B);
    const __nv_bfloat16 *Xg = static_cast<const __nv_bfloat16 *>(a.x);
    const __nv_bfloat16 *Zg = static_cast<const __nv_bfloat16 *>(a.z);
    __nv_bfloat16 *Og = static_cast<__nv_bfloat16 *>(a.out);
    double *lam = reinterpret_cast<double *>(sm + kOffLam);   // first double, then (hi, lo)
    float2 *lam2 = reinterpret_cast<float2 *>(sm + kOffLam);
    float *sdt = reinterpret_cast<float *>(sm + kOffDt);
    float *spt = reinterpret_cast<float *>(sm + kOffPt);
    float *swl = reinterpret_cast<float *>(sm + kOffWl);
    double *stot = reinterpret_cast<double *>(sm + kOffTot);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kOffBar);
    uint32_t *tptr = reinterpret_cast<uint32_t *>(sm + kOffTptr);

    if (warp == 0)
        tmem_alloc(tptr, kCols);
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tptr;
    const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16);   // this warp's lanes

    // ---- the chunk's C and B rows, then its x rows, into shared memory (two commit
    // groups, waited for together); rows past the chunk are zero
    const int nchunks = (L + kL - 1) / kL;
    const int xch = rows / 8;                 // 16-byte chunks of a token's x row
    auto load_cb = [&](int c) {
        const int t0 = c * kL, nt = min(kL, L - t0);
        for (int k = tid; k < kL * 16; k += kThr) {
            const int t = k >> 4, ch = k & 15;
            uint8_t *dc = sm + kOffC + sw128_off(t, ch, kBlkM);
            uint8_t *db = sm + kOffB + sw128_off(t, ch, kBlkM);
            if (t < nt) {
                const int64_t off = (((int64_t)b * T + t0 + t) * G + g) * kNS + ch * 8;
                cp_async16(dc, Cg + off);
                cp_async16(db, Bg + off);
            } else {
                zero16(dc);
                zero16(db);
            }
        }
        cp_async_commit();
    };
    auto load_x = [&](int c) {
        const int t0 = c * kL, nt = min(kL, L - t0);
        for (int k = tid; k < kL * 8; k += kThr) {
            const int t = k >> 3, ch = k & 7;
            uint8_t *dx = sm + kOffXL + t * 128 + ch * 16;
            if (t < nt && ch < xch)
                cp_async16(dx, Xg + (((int64_t)b * T + t0 + t) * H + h) * Dm + row0 + ch * 8);
            else
                zero16(dx);
        }
        cp_async_commit();
    };

    // ---- the state: thread (n = r, half) holds s[d][n] for d = 32 half .. + 31
    S *sbase = static_cast<S *>(a.state) + (int64_t)slot * a.slot_stride +
               ((int64_t)h * Dm + row0) * kNS;
    float st[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int d = 32 * half + j;
        st[j] = d < rows ? ld_f32(sbase, StateCode<S>::v, (int64_t)d * kNS + r) : 0.f;
    }
    // its three pieces, the B operand of D1 (rows d, K = n)
    auto put_state = [&]() {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int d = 32 * half + j;
            __nv_bfloat16 p[kPS];
            split1<kPS>(st[j], p);
            uint8_t *dst = sm + kOffS + (r & 7) * 2;
#pragma unroll
            for (int k = 0; k < kPS; ++k)
                *reinterpret_cast<__nv_bfloat16 *>(dst + sw128_off(k * kDT + d, r >> 3, kPS * kBlkN)) =
                    p[k];
        }
    };
    put_state();
    load_cb(0);
    load_x(0);

    constexpr uint32_t kI64 = idesc_bf16_f32(kL, 64);
    constexpr uint32_t kI192 = idesc_bf16_f32(kL, 3 * kDT);
    constexpr uint32_t kI128 = idesc_bf16_f32(kL, 128);
    const uint32_t base = smem_u32(sm);
    uint32_t ph0 = 0, ph1 = 0;
    int pending = 0;                      // an MMA batch given up on: 1 (D1, D2) or 2 (D3, D4)
    bool complete = true;

    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * kL, nt = min(kL, L - t0);
        // ---- token scalars: dt_eff, the stash's dA and dt, Lambda (prefix sums, double)
        if (tid < kL) {
            float dte = 0.f;
            double l = 0.0;
            if (tid < nt) {
                const int64_t bth = ((int64_t)b * T + t0 + tid) * H + h;
                dte = effective_dt(a.dt[bth], a.dt_bias, h, a.softplus);
                if (write_head) {
                    pa.st_dA[bth] = expf(Ah * dte);
                    pa.st_dt[bth] = dte;
                }
                l = (double)Ah * (double)dte * kLog2e;
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double v = __shfl_up_sync(0xffffffffu, l, o);
                if (lane >= o)
                    l += v;
            }
            sdt[tid] = dte;
            lam[tid] = l;                     // within the warp; warp offsets added below
            if (lane == 31)
                stot[warp] = l;
        }
        cp_async_wait_all();                  // this chunk's C, B and x rows
        fence_async_smem();                   // ... and the state pieces, for the MMAs
        __syncthreads();
        double lfull = 0.0;
        if (tid < kL) {
            double off = 0.0;
            for (int w = 0; w < warp; ++w)
                off += stot[w];
            lfull = lam[tid] + off;
        }
        __syncthreads();                      // every warp total read
        if (tid < kL) {                       // Lambda_t as hi + lo, hi = fp32(Lambda_t)
            const float hi = (float)lfull;
            lam2[tid] = make_float2(hi, (float)(lfull - (double)hi));
        }
        __syncthreads();                      // Lambda complete

        // ---- phase 1: D1 = C s^T, D2 = C B^T (one thread), while the others copy the x
        // rows out of their landing buffer and build B^T, X^T, the per-token factors and
        // the stash's B
        if (tid == 0 && !fault_tx(kFaultPrefill, -1, c)) {
            tc_fence_after();
            uint32_t acc = 0;
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)                   // the pieces stacked
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    tc_mma_bf16(tmem + kD1, desc_k_sw128(base + kOffC + kb * kBlkM + kk * 32),
                                desc_k_sw128(base + kOffS + kb * (kPS * kBlkN) + kk * 32), kI192,
                                acc);
                    acc = 1;
                }
            acc = 0;
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    tc_mma_bf16(tmem + kD2, desc_k_sw128(base + kOffC + kb * kBlkM + kk * 32),
                                desc_k_sw128(base + kOffB + kb * kBlkM + kk * 32), kI128, acc);
                    acc = 1;
                }
            tc_commit(bar);
        }
        {   // the x rows from their landing buffer to the epilogue's buffer, the 16-byte
            // chunks of row t XOR-swizzled by t % 8: the epilogue's lanes read the same
            // chunk of consecutive rows, which then fall on different bank groups
            const uint4 *src = reinterpret_cast<const uint4 *>(sm + kOffXL);
            uint4 *dst = reinterpret_cast<uint4 *>(sm + kOffX);
#pragma unroll
            for (int k = 0; k < kL * 8 / kThr; ++k) {
                const int e = tid + kThr * k, t = e >> 3;
                dst[t * 8 + ((e & 7) ^ (t & 7))] = src[e];
            }
        }
        {   // B^T: one 8 x 8 block per thread. Within each group of 8 lanes the blocks run
            // along a diagonal (n-blocks a, m-blocks a + s), so that both the reads (rows
            // 8 mb + i, chunk nb) and the writes (rows 8 nb + j, chunk mb) of the 8 lanes
            // fall on 8 different 16-byte bank groups of the swizzled layouts
            const int a8 = tid & 7, s8 = (tid >> 3) & 7, mh = (tid >> 6) & 1, nh = tid >> 7;
            const int nb = 8 * nh + a8, mb = 8 * mh + ((a8 + s8) & 7);
            uint4 in[8], out[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                in[i] = *reinterpret_cast<const uint4 *>(sm + kOffB + sw128_off(8 * mb + i, nb, kBlkM));
            transpose8(in, out);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(sm + kOffBT + sw128_off(8 * nb + j, mb, kBlkM)) = out[j];
        }
        if (tid < 128) {   // X^T: 16 token blocks x 8 dim blocks, on diagonals as above
            const int db = tid & 7, tb = 8 * (tid >> 6) + ((db + (tid >> 3)) & 7);
            uint4 in[8], out[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                in[i] = *reinterpret_cast<const uint4 *>(sm + kOffXL + (8 * tb + i) * 128 +
                                                         db * 16);
            transpose8(in, out);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(sm + kOffXT + sw128_off(8 * db + j, tb, kBlkN)) = out[j];
        } else {           // e^{Lambda_t} and w(last, m) dt_m of every token
            const int t = tid - 128;
            const float2 lt = lam2[t], ll = lam2[nt - 1];
            spt[t] = t < nt ? pow2(lt.x + lt.y) : 0.f;
            swl[t] = t < nt ? pow2((ll.x - lt.x) + (ll.y - lt.y)) * sdt[t] : 0.f;
        }
        if (write_group) {   // the stash's B: the chunk's B rows widened
            for (int k = tid; k < nt * 16; k += kThr) {
                const int m = k >> 4, ch = k & 15;
                float f[8];
                Vec16<__nv_bfloat16>::unpack(
                    *reinterpret_cast<const uint4 *>(sm + kOffB + sw128_off(m, ch, kBlkM)), f);
                float *dst = pa.st_B + (((int64_t)b * T + t0 + m) * G + g) * kNS + ch * 8;
                *reinterpret_cast<float4 *>(dst) = make_float4(f[0], f[1], f[2], f[3]);
                *reinterpret_cast<float4 *>(dst + 4) = make_float4(f[4], f[5], f[6], f[7]);
            }
        }
        {
            const bool ok = mbar_wait(bar, ph0);
            if (__syncthreads_or(!ok)) {      // D1 and D2 never completed: give up
                if (tid == 0 && a.err)
                    atomicOr(a.err, SSU_FLAG_TIMEOUT);
                pending = 1;
                complete = false;
                break;
            }
            ph0 ^= 1u;
        }
        tc_fence_after();

        // ---- phase 2: G from D2 (over C and B) and (w dt X)^T (over the state pieces)
        {   // thread (t = r, half): columns m = 64 half .. + 63 of row t. A warp whose 32
            // rows all lie above those columns (or past the chunk) only writes zeros.
            const int t = r;
            const bool zero = 32 * quarter + 31 < 64 * half || 32 * quarter >= nt;
            if (zero) {
#pragma unroll
                for (int jc = 0; jc < 8; ++jc) {
                    const int o = sw128_off(t, 8 * half + jc, kBlkM);
#pragma unroll
                    for (int k = 0; k < kPG; ++k)
                        zero16(sm + kOffG + k * kPieceG + o);
                }
            } else {
                float cbv[2][32];
                tmem_ld32(tl + kD2 + 64 * half, cbv[0]);
                tmem_ld32(tl + kD2 + 64 * half + 32, cbv[1]);
                const float2 lt = lam2[t];
#pragma unroll
                for (int jc = 0; jc < 8; ++jc) {
                    float gv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int m = 64 * half + 8 * jc + e;
                        const float2 lm = lam2[m];
                        gv[e] = (m <= t && t < nt)
                                    ? cbv[jc >> 2][8 * (jc & 3) + e] *
                                          (pow2((lt.x - lm.x) + (lt.y - lm.y)) * sdt[m])
                                    : 0.f;
                    }
                    uint4 p[kPG];
                    split8<kPG>(gv, p);
                    const int o = sw128_off(t, 8 * half + jc, kBlkM);
#pragma unroll
                    for (int k = 0; k < kPG; ++k)
                        *reinterpret_cast<uint4 *>(sm + kOffG + k * kPieceG + o) = p[k];
                }
            }
        }
        for (int k = tid; k < kDT * 16; k += kThr) {   // (d, 8 tokens) per task
            const int d = k >> 4, ch = k & 15;
            const int o = sw128_off(d, ch, kBlkN);
            float xv[8], v[8];
            Vec16<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4 *>(sm + kOffXT + o), xv);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                v[e] = swl[8 * ch + e] * xv[e];
            uint4 p[kPW];
            split8<kPW>(v, p);
#pragma unroll
            for (int q = 0; q < kPW; ++q)
                *reinterpret_cast<uint4 *>(sm + kOffW + sw128_off(q * kDT + d, ch, kPW * kBlkN)) = p[q];
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- phase 3: D3 = G X, D4 = B^T (w dt X) (one thread)
        if (tid == 0) {
            tc_fence_after();
            uint32_t acc = 0;
#pragma unroll
            for (int p = kPG - 1; p >= 0; --p)
#pragma unroll
                for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        tc_mma_bf16(tmem + kD3,
                                    desc_k_sw128(base + kOffG + p * kPieceG + kb * kBlkM + kk * 32),
                                    desc_k_sw128(base + kOffXT + kb * kBlkN + kk * 32), kI64, acc);
                        acc = 1;
                    }
            acc = 0;
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)                   // the pieces stacked
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    tc_mma_bf16(tmem + kD4, desc_k_sw128(base + kOffBT + kb * kBlkM + kk * 32),
                                desc_k_sw128(base + kOffW + kb * (kPW * kBlkN) + kk * 32), kI192,
                                acc);
                    acc = 1;
                }
            tc_commit(bar + 1);
        }
        // this thread's z values (token r, dims 32 half .. + 31) while the products run
        uint4 zr[4];
        {
            const int64_t xi = (((int64_t)b * T + t0 + r) * H + h) * Dm + row0 + 32 * half;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                zr[q] = (Zg && r < nt && 32 * half + 8 * q < rows)
                            ? *reinterpret_cast<const uint4 *>(Zg + xi + 8 * q)
                            : make_uint4(0u, 0u, 0u, 0u);
        }
        {
            const bool ok = mbar_wait(bar + 1, ph1);
            if (__syncthreads_or(!ok)) {      // D3 and D4 never completed: give up
                if (tid == 0 && a.err)
                    atomicOr(a.err, SSU_FLAG_TIMEOUT);
                pending = 2;
                complete = false;
                break;
            }
            ph1 ^= 1u;
        }
        tc_fence_after();
        if (c + 1 < nchunks) {                // C, B and G (the x landing buffer) are free
            load_cb(c + 1);
            load_x(c + 1);
        }

        // ---- phase 4: outputs of token t = r, dims 32 half .. + 31
        {
            float d1[32], d3[32];
            tmem_ld32(tl + kD1 + 2 * kDT + 32 * half, d1);          // pieces, smallest first
#pragma unroll
            for (int p = kPS - 2; p >= 0; --p) {
                float dp[32];
                tmem_ld32(tl + kD1 + p * kDT + 32 * half, dp);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    d1[j] += dp[j];
            }
            tmem_ld32(tl + kD3 + 32 * half, d3);
            const int t = r;
            if (t < nt) {
                const int64_t xi = (((int64_t)b * T + t0 + t) * H + h) * Dm + row0 + 32 * half;
                const float pt = spt[t];
                float xv[32], y[32];
                const uint8_t *xrow = sm + kOffX + t * 128;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    Vec16<__nv_bfloat16>::unpack(
                        *reinterpret_cast<const uint4 *>(xrow + (((4 * half + q) ^ (t & 7)) << 4)),
                        xv + 8 * q);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    y[j] = fmaf(pt, d1[j], d3[j]) + Dh * xv[j];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (32 * half + 8 * q >= rows)
                        break;
                    if (Zg) {
                        float zf[8];
                        Vec16<__nv_bfloat16>::unpack(zr[q], zf);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            y[8 * q + e] *= __fdividef(zf[e], 1.f + __expf(-zf[e]));
                    }
                    float yy[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        yy[e] = y[8 * q + e];
                    *reinterpret_cast<uint4 *>(Og + xi + 8 * q) = Vec16<__nv_bfloat16>::pack(yy);
                    if (stash) {
                        float *u = pa.st_U + xi + 8 * q;
                        *reinterpret_cast<float4 *>(u) =
                            make_float4(xv[8 * q], xv[8 * q + 1], xv[8 * q + 2], xv[8 * q + 3]);
                        *reinterpret_cast<float4 *>(u + 4) =
                            make_float4(xv[8 * q + 4], xv[8 * q + 5], xv[8 * q + 6], xv[8 * q + 7]);
                    }
                }
            }
        }
        // ---- the state: s[d][n] = e^{Lambda_last} s[d][n] + D4[n][d], then its pieces
        {
            float d4[32];
            tmem_ld32(tl + kD4 + 2 * kDT + 32 * half, d4);          // pieces, smallest first
#pragma unroll
            for (int p = kPW - 2; p >= 0; --p) {
                float dp[32];
                tmem_ld32(tl + kD4 + p * kDT + 32 * half, dp);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    d4[j] += dp[j];
            }
            const float pl = spt[nt - 1];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                st[j] = fmaf(pl, st[j], d4[j]);
            if (c + 1 < nchunks)
                put_state();
        }
        tc_fence_before();
        fence_async_smem();
        __syncthreads();                      // this chunk's x rows and accumulators are read
    }

    // ---- the final state, once (the stash mode leaves the committed state read-only)
    if (complete && !stash) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int d = 32 * half + j;
            if (d < rows)
                st_f32(sbase, StateCode<S>::v, (int64_t)d * kNS + r, st[j]);
        }
    }
    // After a give-up, the MMA batch it gave up on is waited for once more (bounded)
    // before the tensor memory is released; should that wait run out too (never
    // expected), those MMAs may still write the released columns.
    if (pending == 1)
        mbar_wait(bar, ph0);
    else if (pending == 2)
        mbar_wait(bar + 1, ph1);
    cp_async_wait_all();                      // no copy outlives the CTA
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        tmem_dealloc(tmem, kCols);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

template <typename S>
int launch_s(const PrefillArgs &a, cudaStream_t stream)
{
    const int dtiles = (a.d.Dm + kDT - 1) / kDT;
    const int64_t grid = (int64_t)a.d.active * a.d.H * dtiles;
    if (grid == 0 || a.T == 0)
        return SSU_OK;
    if (grid > 0x7fffffffLL)
        return SSU_ERR_SHAPE;
    const KernelFacts *f = kernel_facts<ssu_prefill_tc_kernel<S>>(kThr, kSmem);
    if (!f || f->status != SSU_OK)
        return SSU_ERR_CUDA;
    return launch_kernel(ssu_prefill_tc_kernel<S>, (unsigned)grid, kThr, kSmem, stream, a,
                         dtiles);
}

}  // namespace

#ifdef SSU_WAIT_TEST
SSU_WAIT_FAULT_SETTER(wait_fault_set_prefill_tc)
#endif

// The chunked tensor-core form when it applies (bf16 x, z, B and C; dstate 128; dim a
// multiple of 8; 16-byte aligned rows of x, z, out and the stash's U); -1 otherwise.
int launch_prefill_tc(const PrefillArgs &a, int state_dtype, cudaStream_t s)
{
    const DecodeArgs &d = a.d;
    if (d.N != kNS || d.x_dtype != SSU_BF16 || d.bc_dtype != SSU_BF16 || d.Dm % 8 != 0)
        return -1;
    if (!aligned16(d.x) || !aligned16(d.out) || !aligned16(d.B) || !aligned16(d.C) ||
        (d.z && !aligned16(d.z)) || (a.st_U && !aligned16(a.st_U)) ||
        (a.st_B && !aligned16(a.st_B)))
        return -1;
    switch (state_dtype) {
    case SSU_F32: return launch_s<float>(a, s);
    case SSU_F16: return launch_s<__half>(a, s);
    case SSU_BF16: return launch_s<__nv_bfloat16>(a, s);
    default: return SSU_ERR_DTYPE;
    }
}

}  // namespace ssu
