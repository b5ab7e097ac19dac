// ssu_ddtree.cu -- tree verify: the output of every node of a draft tree, each from the
// committed state along its own ancestor path, in one launch.
//
// Selective State Update page (TensorRT-Edge-LLM C++ API),
// mamba_ssm::invokeSelectiveStateUpdateDDTree: the committed state stays read-only; for
// every verify node the recurrence runs from the committed state over the node's
// ancestor path in root-to-node order, the node's output is taken there, and the node's
// own (dA, x, B, dt) tuple goes to the replay stash for the accepted-path commit. Trees
// hold at most 128 nodes.
//
// Walking every path separately would cost one full state update per path node. The
// kernel unrolls the recurrence along the path j_0 .. j_k = i instead:
//     s_i = W_i * s0 + sum_m w_im * dt_jm * x_jm * B_jm,
//     w_im = product of dA_jl over l > m,   W_i = product of dA over the whole path,
// so that with a_i = s0 . C_i (one dot product over dstate per dim row)
//     out_i = W_i * a_i + sum_m w_im * dt_jm * (C_i . B_jm) * x_jm + D * x_i.
// The only dense work is a_i, dim x dstate multiply-adds per node and head (one decode
// step without its state write); the path sums cost (path length) x (dim + dstate). No
// node's state is ever formed and nothing is written to the pool.
//
// Work items are (row, head, 64-row dim tile), row-major. A persistent CTA of 8 warps
// takes a contiguous range of items, so consecutive items share their row's tree and its
// C . B products, built once per (row, group) in shared memory:
//   * parents of the row, each node's path checked (exactly depth parent steps, then
//     parent -1; otherwise the node is malformed: outputs 0, SSU_FLAG_TREE);
//   * C of every node widened to fp32 (rows padded against bank conflicts);
//   * for every node i and every node j_m on its path: j_m and cb = C_i . B_jm.
// Per item, the path coefficients w_im * dt_jm * cb and W_i are formed once per node;
// a lane holds two dim rows of the committed state over one column group (64 columns at
// dstate 128) in registers and accumulates a_i with packed FP32 FMAs against broadcast
// shared loads of C_i; the column groups' partial sums meet in shared memory, and the
// epilogue adds the path sums and writes the outputs.
#include "ssu_common.cuh"

namespace ssu {
namespace {

constexpr int kThreads = 256;      // 8 warps, one CTA per SM
constexpr int kTile = 64;          // dim rows per work item, two per lane
constexpr int kMaxNodes = 128;     // the verify budget
constexpr int kChunk = 16;         // nodes whose a_i are formed between two barriers

template <int N> struct TGeo {
    static constexpr int CH = N > 64 ? N / 64 : 1;    // column groups
    static constexpr int K = N / CH;                  // state columns per lane
    static constexpr int NG = (kThreads / 32) / CH;   // node groups
    static constexpr int NPG = kChunk / NG;           // nodes per group and chunk
    static constexpr int CP = N + 4;                  // padded fp32 row of C (floats)
    static_assert(K % 4 == 0 && NPG >= 1 && NG * NPG == kChunk, "tree geometry");
};

// Shared-memory layout (byte offsets, 16-byte aligned). E = T (T + 1) / 2 bounds the
// number of (node, path node) pairs.
struct TLayout {
    int cf, xs, cb, coef, pj, part, par, cnt, off, da, dtv, wt, total;
    __host__ __device__ static int up16(int v) { return (v + 15) & ~15; }
    __host__ __device__ TLayout(int T, int N, int ch, int es_x)
    {
        const int E = T * (T + 1) / 2;
        cf = 0;
        xs = cf + up16(T * (N + 4) * 4);
        cb = xs + up16(T * kTile * es_x);
        coef = cb + up16(E * 4);
        pj = coef + up16(E * 4);
        part = pj + up16(E * 2);
        par = part + ch * kChunk * kTile * 4;
        cnt = par + up16(T * 4);
        off = cnt + up16(T * 4);
        da = off + up16(T * 4);
        dtv = da + up16(T * 4);
        wt = dtv + up16(T * 4);
        total = wt + up16(T * 4);
    }
};

// C_i . B_j over dstate: C_i from shared memory (fp32), B_j from global memory (16-byte
// rows of the input type).
template <int N>
__device__ __forceinline__ float dot_cb(const float *ci, const void *B, int dtype,
                                        int64_t base)
{
    float s0 = 0.f, s1 = 0.f;
    if (dtype == SSU_F32) {
        const float4 *bp = reinterpret_cast<const float4 *>(static_cast<const float *>(B) + base);
#pragma unroll 4
        for (int q = 0; q < N / 4; ++q) {
            const float4 bv = __ldg(bp + q);
            const float4 cv = *reinterpret_cast<const float4 *>(ci + 4 * q);
            s0 = fmaf(cv.x, bv.x, s0);
            s1 = fmaf(cv.y, bv.y, s1);
            s0 = fmaf(cv.z, bv.z, s0);
            s1 = fmaf(cv.w, bv.w, s1);
        }
    } else {
        const uint4 *bp =
            reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(B) + base);
#pragma unroll 2
        for (int q = 0; q < N / 8; ++q) {
            const uint4 raw = __ldg(bp + q);
            float f[8];
            if (dtype == SSU_BF16)
                Vec16<__nv_bfloat16>::unpack(raw, f);
            else
                Vec16<__half>::unpack(raw, f);
            const float4 c0 = *reinterpret_cast<const float4 *>(ci + 8 * q);
            const float4 c1 = *reinterpret_cast<const float4 *>(ci + 8 * q + 4);
            s0 = fmaf(c0.x, f[0], s0);
            s1 = fmaf(c0.y, f[1], s1);
            s0 = fmaf(c0.z, f[2], s0);
            s1 = fmaf(c0.w, f[3], s1);
            s0 = fmaf(c1.x, f[4], s0);
            s1 = fmaf(c1.y, f[5], s1);
            s0 = fmaf(c1.z, f[6], s0);
            s1 = fmaf(c1.w, f[7], s1);
        }
    }
    return s0 + s1;
}

// Element e of the x tile held in shared memory in its input type.
__device__ __forceinline__ float xs_at(const uint8_t *xs, int x_dtype, int e)
{
    if (x_dtype == SSU_F32)
        return reinterpret_cast<const float *>(xs)[e];
    return bits_f32(reinterpret_cast<const uint16_t *>(xs)[e], x_dtype);
}

// Shared state of one (row, group): parents, path checks, C, path nodes and C . B.
template <int N>
__device__ void stage_row(const TreeArgs &ta, const TLayout &lay, uint8_t *sm, int b, int g,
                          bool reporter)
{
    using Gm = TGeo<N>;
    const DecodeArgs &a = ta.d;
    const int T = ta.T, G = a.G, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *Cf = reinterpret_cast<float *>(sm + lay.cf);
    float *cb = reinterpret_cast<float *>(sm + lay.cb);
    uint16_t *pj = reinterpret_cast<uint16_t *>(sm + lay.pj);
    int *par = reinterpret_cast<int *>(sm + lay.par);
    int *cnt = reinterpret_cast<int *>(sm + lay.cnt);
    int *off = reinterpret_cast<int *>(sm + lay.off);

    for (int i = tid; i < T; i += kThreads)
        par[i] = ta.parents[(int64_t)b * T + i];
    for (int e = tid; e < T * N; e += kThreads) {
        const int i = e / N, n = e % N;
        Cf[i * Gm::CP + n] = ld_f32(a.C, a.bc_dtype, (((int64_t)b * T + i) * G + g) * N + n);
    }
    __syncthreads();
    // every node's walk: exactly depth parent steps inside [0, T), then parent -1
    for (int i = tid; i < T; i += kThreads) {
        const int depth = ta.depths[(int64_t)b * T + i];
        bool ok = depth >= 0 && depth < kMaxNodes;
        int j = i;
        for (int k = 0; ok && k < depth; ++k) {
            j = par[j];
            ok = j >= 0 && j < T;
        }
        ok = ok && par[j] == -1;
        cnt[i] = ok ? depth + 1 : 0;
        if (!ok && reporter && a.err)
            atomicOr(a.err, SSU_FLAG_TREE);
    }
    __syncthreads();
    if (warp == 0) {                     // exclusive prefix sum of the path lengths
        int carry = 0;
        for (int base = 0; base < T; base += 32) {
            const int i = base + lane;
            const int v = i < T ? cnt[i] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += t;
            }
            if (i < T)
                off[i] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    __syncthreads();
    // path nodes and C_i . B_j: two threads per node, alternate path entries
    for (int t = tid; t < 2 * T; t += kThreads) {
        const int i = t >> 1, p = t & 1, c = cnt[i], o = off[i];
        int j = i;
        for (int k = 0; k < c; ++k) {
            if ((k & 1) == p) {
                pj[o + k] = static_cast<uint16_t>(j);
                cb[o + k] = dot_cb<N>(Cf + i * Gm::CP, a.B, a.bc_dtype,
                                      (((int64_t)b * T + j) * G + g) * N);
            }
            j = par[j];
        }
    }
}

// Per-item values: dt_eff and dA of every node for head h (and their stash entries), the
// x tile (and the U stash), the B stash once per (row, group).
__device__ void stage_item(const TreeArgs &ta, const TLayout &lay, uint8_t *sm, int b, int h,
                           int g, int row0, int rows, int dtile)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, G = a.G, Dm = a.Dm, N = a.N, tid = threadIdx.x;
    const int es_x = a.x_dtype == SSU_F32 ? 4 : 2;
    uint8_t *Xs = sm + lay.xs;
    float *sdA = reinterpret_cast<float *>(sm + lay.da);
    float *sdt = reinterpret_cast<float *>(sm + lay.dtv);
    const float Ah = a.A[h];
    for (int i = tid; i < T; i += kThreads) {
        const int64_t bi = (int64_t)b * T + i;
        const float dte = effective_dt(a.dt[bi * H + h], a.dt_bias, h, a.softplus);
        const float dA = expf(Ah * dte);
        sdA[i] = dA;
        sdt[i] = dte;
        if (dtile == 0) {
            ta.st_dA[bi * H + h] = dA;
            ta.st_dt[bi * H + h] = dte;
        }
    }
    for (int e = tid; e < T * kTile; e += kThreads) {
        const int i = e / kTile, d = e % kTile;
        uint32_t v = 0;
        if (d < rows) {
            const int64_t xi = (((int64_t)b * T + i) * H + h) * Dm + row0 + d;
            v = ld_bits(a.x, a.x_dtype, xi);
            ta.st_U[xi] = bits_f32(v, a.x_dtype);
        }
        if (es_x == 4)
            reinterpret_cast<uint32_t *>(Xs)[e] = v;
        else
            reinterpret_cast<uint16_t *>(Xs)[e] = static_cast<uint16_t>(v);
    }
    if (dtile == 0 && h % (H / G) == 0) {
        for (int e = tid; e < T * N; e += kThreads) {
            const int64_t bi = ((int64_t)b * T + e / N) * G + g;
            ta.st_B[bi * N + e % N] = ld_f32(a.B, a.bc_dtype, bi * N + e % N);
        }
    }
}

// Path coefficients of head h: coef[o_i + m] = w_im * dt_jm * cb[o_i + m], W_i.
__device__ void path_coefs(const TLayout &lay, uint8_t *sm, int T)
{
    const float *cb = reinterpret_cast<const float *>(sm + lay.cb);
    float *coef = reinterpret_cast<float *>(sm + lay.coef);
    const uint16_t *pj = reinterpret_cast<const uint16_t *>(sm + lay.pj);
    const int *cnt = reinterpret_cast<const int *>(sm + lay.cnt);
    const int *off = reinterpret_cast<const int *>(sm + lay.off);
    const float *sdA = reinterpret_cast<const float *>(sm + lay.da);
    const float *sdt = reinterpret_cast<const float *>(sm + lay.dtv);
    float *wt = reinterpret_cast<float *>(sm + lay.wt);
    for (int i = threadIdx.x; i < T; i += kThreads) {
        const int c = cnt[i], o = off[i];
        float w = 1.f;
        for (int k = 0; k < c; ++k) {
            const int j = pj[o + k];
            coef[o + k] = w * sdt[j] * cb[o + k];
            w *= sdA[j];
        }
        wt[i] = w;
    }
}

template <typename S, int N>
__global__ void __launch_bounds__(kThreads, 1)
ssu_ddtree_kernel(const __grid_constant__ TreeArgs ta, const int dtiles, const int64_t nitems)
{
    using Gm = TGeo<N>;
    extern __shared__ __align__(16) uint8_t sm[];
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, Dm = a.Dm, hpg = H / a.G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ch = warp % Gm::CH, ng = warp / Gm::CH;
    const int es_x = a.x_dtype == SSU_F32 ? 4 : 2;
    const TLayout lay(T, N, Gm::CH, es_x);
    const float *Cf = reinterpret_cast<const float *>(sm + lay.cf);
    const uint8_t *Xs = sm + lay.xs;
    const float *coef = reinterpret_cast<const float *>(sm + lay.coef);
    const uint16_t *pj = reinterpret_cast<const uint16_t *>(sm + lay.pj);
    float *part = reinterpret_cast<float *>(sm + lay.part);
    const int *cnt = reinterpret_cast<const int *>(sm + lay.cnt);
    const int *off = reinterpret_cast<const int *>(sm + lay.off);
    const float *wt = reinterpret_cast<const float *>(sm + lay.wt);

    const int64_t first = nitems * blockIdx.x / gridDim.x;
    const int64_t last = nitems * (blockIdx.x + 1) / gridDim.x;
    int cur_b = -1, cur_g = -1;
    for (int64_t it = first; it < last; ++it) {
        const int dtile = (int)(it % dtiles);
        const int h = (int)((it / dtiles) % H);
        const int b = (int)(it / ((int64_t)dtiles * H));
        const int g = h / hpg;
        const int row0 = dtile * kTile;
        const int rows = min(kTile, Dm - row0);
        const bool reporter = h == 0 && dtile == 0;
        const int slot = a.idx ? a.idx[b] : b;
        if (slot < 0) {                  // padding row: zero outputs at every node
            for (int e = tid; e < T * rows; e += kThreads) {
                const int i = e / rows, d = e % rows;
                st_f32(a.out, a.x_dtype, (((int64_t)b * T + i) * H + h) * Dm + row0 + d, 0.f);
            }
            continue;
        }
        if (slot >= a.P) {
            if (reporter && tid == 0 && a.err)
                atomicOr(a.err, SSU_FLAG_INDEX_RANGE);
            continue;
        }
        __syncthreads();                 // shared memory of the previous item is free
        if (b != cur_b || g != cur_g) {
            stage_row<N>(ta, lay, sm, b, g, reporter);
            cur_b = b;
            cur_g = g;
        }
        stage_item(ta, lay, sm, b, h, g, row0, rows, dtile);

        // the lane's two dim rows of the committed state, one column group
        const S *base = static_cast<const S *>(a.state) + (int64_t)slot * a.slot_stride +
                        (int64_t)h * Dm * N + ch * Gm::K;
        float2 s[2][Gm::K / 2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int d = lane + 32 * r;
#pragma unroll
            for (int q = 0; q < Gm::K / 4; ++q) {
                const float4 v = d < rows ? Quad<S>::load(base + (int64_t)(row0 + d) * N + 4 * q)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                s[r][2 * q] = make_float2(v.x, v.y);
                s[r][2 * q + 1] = make_float2(v.z, v.w);
            }
        }
        __syncthreads();                 // sdA, sdt, x tile (and the row's tables) ready
        path_coefs(lay, sm, T);
        const float Dh = a.D ? a.D[h] : 0.f;

        const int nchunks = (T + kChunk - 1) / kChunk;
        for (int c = 0; c < nchunks; ++c) {
            // ---- a_i over this warp's column group for its NPG nodes of the chunk
            const int n0 = c * kChunk + ng * Gm::NPG;
            const float *crow[Gm::NPG];
#pragma unroll
            for (int nd = 0; nd < Gm::NPG; ++nd)
                crow[nd] = Cf + (n0 + nd < T ? n0 + nd : 0) * Gm::CP + ch * Gm::K;
            float2 acc[Gm::NPG][2];
#pragma unroll
            for (int nd = 0; nd < Gm::NPG; ++nd)
                acc[nd][0] = acc[nd][1] = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < Gm::K / 4; ++q) {
#pragma unroll
                for (int nd = 0; nd < Gm::NPG; ++nd) {
                    const float4 cv = *reinterpret_cast<const float4 *>(crow[nd] + 4 * q);
                    const float2 lo = make_float2(cv.x, cv.y), hi = make_float2(cv.z, cv.w);
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        acc[nd][r] = __ffma2_rn(s[r][2 * q], lo, acc[nd][r]);
                        acc[nd][r] = __ffma2_rn(s[r][2 * q + 1], hi, acc[nd][r]);
                    }
                }
            }
#pragma unroll
            for (int nd = 0; nd < Gm::NPG; ++nd)
#pragma unroll
                for (int r = 0; r < 2; ++r)
                    part[(ch * kChunk + ng * Gm::NPG + nd) * kTile + lane + 32 * r] =
                        acc[nd][r].x + acc[nd][r].y;
            __syncthreads();                 // partial sums (and path coefficients) ready

            // ---- epilogue: out_i = W_i a_i + sum over the path + D x_i
            for (int e = tid; e < kChunk * kTile; e += kThreads) {
                const int n = e / kTile, d = e % kTile, i = c * kChunk + n;
                if (i >= T || d >= rows)
                    continue;
                float av = 0.f;
#pragma unroll
                for (int q = 0; q < Gm::CH; ++q)
                    av += part[(q * kChunk + n) * kTile + d];
                float y = 0.f;
                const int cn = cnt[i];
                if (cn > 0) {
                    const int o = off[i];
                    float p0 = 0.f, p1 = 0.f;
                    int k = 0;
                    for (; k + 1 < cn; k += 2) {
                        p0 = fmaf(coef[o + k], xs_at(Xs, a.x_dtype, pj[o + k] * kTile + d), p0);
                        p1 = fmaf(coef[o + k + 1],
                                  xs_at(Xs, a.x_dtype, pj[o + k + 1] * kTile + d), p1);
                    }
                    if (k < cn)
                        p0 = fmaf(coef[o + k], xs_at(Xs, a.x_dtype, pj[o + k] * kTile + d), p0);
                    y = fmaf(wt[i], av, p0 + p1) + Dh * xs_at(Xs, a.x_dtype, i * kTile + d);
                }
                st_f32(a.out, a.x_dtype, (((int64_t)b * T + i) * H + h) * Dm + row0 + d, y);
            }
            __syncthreads();                 // part is free for the next chunk
        }
    }
}

template <typename S, int N>
int launch_n(const TreeArgs &a, cudaStream_t stream)
{
    using Gm = TGeo<N>;
    const int dtiles = (a.d.Dm + kTile - 1) / kTile;
    const int64_t nitems = (int64_t)a.d.active * a.d.H * dtiles;
    if (nitems == 0 || a.T == 0)
        return SSU_OK;
    const int es_x = a.d.x_dtype == SSU_F32 ? 4 : 2;
    const TLayout lay(a.T, N, Gm::CH, es_x);
    if (lay.total > 227 * 1024)
        return SSU_ERR_UNSUPPORTED;
    static int configured[64], sms[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        dev = 0;
    if (configured[dev] < lay.total) {
        if (cudaFuncSetAttribute(ssu_ddtree_kernel<S, N>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 227 * 1024) != cudaSuccess)
            return SSU_ERR_CUDA;
        configured[dev] = 227 * 1024;
    }
    if (sms[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        sms[dev] = n > 0 ? n : 148;
    }
    const int64_t grid = nitems < sms[dev] ? nitems : sms[dev];
    ssu_ddtree_kernel<S, N><<<(unsigned)grid, kThreads, lay.total, stream>>>(a, dtiles, nitems);
    return SSU_OK;
}

template <typename S>
int launch_s(const TreeArgs &a, cudaStream_t s)
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

int launch_ddtree(const TreeArgs &a, int state_dtype, cudaStream_t s)
{
    switch (state_dtype) {
    case SSU_F32: return launch_s<float>(a, s);
    case SSU_F16: return launch_s<__half>(a, s);
    case SSU_BF16: return launch_s<__nv_bfloat16>(a, s);
    default: return SSU_ERR_DTYPE;
    }
}

}  // namespace ssu
